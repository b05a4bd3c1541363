"""Seeded synthetic video-token workloads for block-sparse Top-p attention.

This module only draws random tensors; it holds none of the method's arithmetic
(no pooling, scoring, softmax, selection or attention). Both the CPU oracle and
the CUDA path consume the tensors it returns.

Structure of the inputs (per the workloads the pages describe: video DiT layers whose
latent frames are rasters of tokens, FVAttn page "AI视频生成的阿喀琉斯之踵" section):

    Q[b,h,t,:] = tau_h * (N_Q + alpha_h * c[frame(t), region(t)])
    K[b,h,t,:] =          N_K + alpha_h * c[frame(t), region(t)]
    V[b,h,t,:] = N_V

with N_* i.i.d. standard normal, frame(t) = t // frame_len, region(t) = (t mod frame_len) //
region_len, and one centroid c ~ N(0, I_d) per (frame, region), shared by Q, K and all heads.
alpha_h and tau_h are per-head draws (or constants). Draw order is fixed: N_Q, N_K, N_V,
centroids, alpha, tau. Generation can run on the CPU or on a CUDA device (torch Philox);
the two give different but individually reproducible values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import torch

__all__ = ["Workload", "WORKLOADS", "get_workload", "make_inputs", "P_SWEEP"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    d: int
    frame_len: int
    region_len: int
    dtype: str                      # "f32" or "bf16"
    alpha: Tuple                    # ("const", a) or ("uniform", lo, hi)
    tau: Optional[Tuple] = None     # None or ("logu", lo, hi)
    seed: int = 0
    p: float = 0.9
    block: int = 64

    @property
    def frames(self) -> int:
        return -(-self.S // self.frame_len)

    @property
    def nb(self) -> int:
        return -(-self.S // self.block)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the layer study. Sizes: tokens per latent frame are given by the
# latent raster (30x52 = 1560, 45x80 = 3600).
WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=2, S=1024, d=64, frame_len=256, region_len=64,
                     dtype="f32", alpha=("const", 2.0), seed=0),
    "single": Workload("single", B=1, H=12, S=8192, d=128, frame_len=1024, region_len=256,
                       dtype="bf16", alpha=("uniform", 0.0, 3.0), seed=1),
    "dit": Workload("dit", B=1, H=40, S=32760, d=128, frame_len=1560, region_len=256,
                    dtype="bf16", alpha=("uniform", 0.0, 3.0), tau=("logu", 0.5, 4.0), seed=2),
    "psweep": Workload("psweep", B=1, H=12, S=32760, d=128, frame_len=1560, region_len=256,
                       dtype="bf16", alpha=("uniform", 0.0, 3.0), seed=3),
    "long": Workload("long", B=1, H=40, S=75600, d=128, frame_len=3600, region_len=256,
                     dtype="bf16", alpha=("uniform", 0.0, 3.0), seed=4),
}

P_SWEEP = (0.5, 0.8, 0.9, 0.95, 0.99, 1.0)


def get_workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.replace(**overrides) if overrides else w


def _torch_dtype(s: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[s]


def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None):
    """Draw (Q, K, V) of shape [B, H, S, d] in w.dtype on `device`, plus the per-head draws.

    Returns a dict with q, k, v (contiguous), alpha [H] and tau [H] (fp32, on the CPU).
    """
    seed = w.seed if seed is None else seed
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    shape = (w.B, w.H, w.S, w.d)
    f32 = torch.float32
    nq = torch.randn(shape, generator=g, device=dev, dtype=f32)
    nk = torch.randn(shape, generator=g, device=dev, dtype=f32)
    v = torch.randn(shape, generator=g, device=dev, dtype=f32)
    regions = -(-w.frame_len // w.region_len)
    cent = torch.randn((w.frames, regions, w.d), generator=g, device=dev, dtype=f32)
    if w.alpha[0] == "const":
        alpha = torch.full((w.H,), float(w.alpha[1]), device=dev, dtype=f32)
    elif w.alpha[0] == "uniform":
        lo, hi = w.alpha[1], w.alpha[2]
        alpha = lo + (hi - lo) * torch.rand((w.H,), generator=g, device=dev, dtype=f32)
    else:
        raise ValueError(w.alpha)
    if w.tau is None:
        tau = torch.ones((w.H,), device=dev, dtype=f32)
    elif w.tau[0] == "logu":
        lo, hi = math.log(w.tau[1]), math.log(w.tau[2])
        tau = torch.exp(lo + (hi - lo) * torch.rand((w.H,), generator=g, device=dev, dtype=f32))
    else:
        raise ValueError(w.tau)

    t = torch.arange(w.S, device=dev)
    fr = t // w.frame_len
    rg = (t % w.frame_len) // w.region_len
    c_tok = cent[fr, rg]                                   # [S, d]
    a = alpha.view(1, w.H, 1, 1)
    struct = a * c_tok.view(1, 1, w.S, w.d)                # [1, H, S, d]
    q = (nq + struct) * tau.view(1, w.H, 1, 1)
    k = nk + struct
    del nq, nk, struct
    dt = _torch_dtype(w.dtype)
    return {
        "q": q.to(dt).contiguous(),
        "k": k.to(dt).contiguous(),
        "v": v.to(dt).contiguous(),
        "alpha": alpha.cpu(),
        "tau": tau.cpu(),
    }
