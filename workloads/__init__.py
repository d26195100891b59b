"""Seeded synthetic inputs for the KDA core.

This module is shared by the CUDA path's tests/bench and by the oracle's tests.
It holds none of the method's arithmetic: it only draws random numbers, in a
fixed order, and rounds them to the input dtype.  Every normalisation,
sigmoid and gate is applied by the library's in-kernel switches on the GPU and,
independently, by the oracle in float64.

Workloads (sizes from the KDA layer geometry Dk = Dv = 128 of Kimi K3):
  tiny_fp32      B=1  H=HV=2   T=64     D=16  C=16  fp32, A_log=0, S0=0, seed 0
  prefill_bf16   B=1  H=HV=16  T=4096   D=128 C=64  bf16, A_log~U(-1,1), S0~N(0,0.02)
  gva_bf16       B=4  H=16 HV=32 T=8192 D=128 C=64  bf16, A_log~U(-1,1), dt_bias~N(0,0.5)
  kcp_bf16       B=1  H=HV=16  T=65536 (8 x 8192) D=128 C=64 bf16, as prefill
  decode_bf16    B=256 H=HV=32 D=128, S~N(0,0.05) fp32, 512 steps, bf16 q/k/v

Draw order: q, k, v, z, beta-logit, A_log, dt_bias, S0 (one torch.Generator per
workload, seeded with the workload index unless stated).  N(0, s) means standard
deviation s.  q, k, v, z and beta-logits are N(0,1) unless a caller overrides
their distribution for an edge case.
"""
from dataclasses import dataclass, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    HV: int
    Dk: int
    Dv: int
    chunk: int
    dtype: str            # "f32" or "bf16": dtype of q, k, v, z, beta and o
    seed: int
    a_log: str = "zero"   # "zero" or "uniform" (U(-1,1) per value head)
    dt_bias_std: Optional[float] = None
    s0_std: Optional[float] = None
    n_seg: int = 1
    steps: int = 0        # decode workloads: consecutive steps

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def token_heads(self) -> int:
        return self.B * self.T * self.HV


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", B=1, T=64, H=2, HV=2, Dk=16, Dv=16, chunk=16,
                          dtype="f32", seed=0),
    "prefill_bf16": Workload("prefill_bf16", B=1, T=4096, H=16, HV=16, Dk=128, Dv=128,
                             chunk=64, dtype="bf16", seed=1, a_log="uniform", s0_std=0.02),
    "gva_bf16": Workload("gva_bf16", B=4, T=8192, H=16, HV=32, Dk=128, Dv=128, chunk=64,
                         dtype="bf16", seed=2, a_log="uniform", dt_bias_std=0.5),
    "kcp_bf16": Workload("kcp_bf16", B=1, T=65536, H=16, HV=16, Dk=128, Dv=128, chunk=64,
                         dtype="bf16", seed=3, a_log="uniform", s0_std=0.02, n_seg=8),
    "decode_bf16": Workload("decode_bf16", B=256, T=1, H=32, HV=32, Dk=128, Dv=128, chunk=1,
                            dtype="bf16", seed=4, s0_std=0.05, steps=512),
}
ORDER = ["tiny_fp32", "prefill_bf16", "gva_bf16", "kcp_bf16", "decode_bf16"]


def workload(name: str, **overrides) -> Workload:
    """A named workload, optionally with fields replaced (e.g. a smaller T)."""
    return replace(WORKLOADS[name], **overrides) if overrides else WORKLOADS[name]


def _normal(gen, shape, std=1.0, mean=0.0, device="cpu"):
    x = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x


def _uniform(gen, shape, lo, hi, device="cpu"):
    x = torch.rand(shape, generator=gen, dtype=torch.float32, device=device)
    return x.mul_(hi - lo).add_(lo)


def chunk_inputs(w: Workload, seed: Optional[int] = None, device="cpu",
                 z_mean: float = 0.0, z_std: float = 1.0):
    """Raw inputs for one chunked forward of workload ``w``.

    Returns a dict of tensors on ``device``:
      q, k [B,T,H,Dk], v [B,T,HV,Dv], g (raw gate input z) [B,T,HV,Dk],
      beta (logit) [B,T,HV]  -- all in w's dtype;
      A_log [HV] fp32, dt_bias [HV,Dk] fp32 or None, S0 [B,HV,Dk,Dv] fp32 or None.
    All three in-kernel switches are meant to be on for these inputs.
    ``z_mean``/``z_std`` shift the gate input (slow- or fast-decay edge cases).
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed if seed is None else seed)
    dt = w.torch_dtype
    B, T, H, HV, Dk, Dv = w.B, w.T, w.H, w.HV, w.Dk, w.Dv
    q = _normal(gen, (B, T, H, Dk), device=device).to(dt)
    k = _normal(gen, (B, T, H, Dk), device=device).to(dt)
    v = _normal(gen, (B, T, HV, Dv), device=device).to(dt)
    z = _normal(gen, (B, T, HV, Dk), std=z_std, mean=z_mean, device=device).to(dt)
    beta = _normal(gen, (B, T, HV), device=device).to(dt)
    if w.a_log == "uniform":
        A_log = _uniform(gen, (HV,), -1.0, 1.0, device=device)
    else:
        A_log = torch.zeros(HV, dtype=torch.float32, device=device)
    dt_bias = (_normal(gen, (HV, Dk), std=w.dt_bias_std, device=device)
               if w.dt_bias_std is not None else None)
    S0 = (_normal(gen, (B, HV, Dk, Dv), std=w.s0_std, device=device)
          if w.s0_std is not None else None)
    return {"q": q, "k": k, "v": v, "g": z, "beta": beta, "A_log": A_log,
            "dt_bias": dt_bias, "S0": S0}


def activated_inputs(w: Workload, seed: Optional[int] = None, device="cpu", g_min=-5.0):
    """Inputs for the switches-off path: values drawn directly in the ranges the
    switches would produce, with no arithmetic of the method applied.

      q, k ~ N(0, 1/Dk) (near-unit norm), v ~ N(0,1),
      g ~ U(g_min, 0) (log-decay), beta ~ U(0,1), S0 as the workload says.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed if seed is None else seed)
    dt = w.torch_dtype
    B, T, H, HV, Dk, Dv = w.B, w.T, w.H, w.HV, w.Dk, w.Dv
    s = 1.0 / (Dk ** 0.5)
    q = _normal(gen, (B, T, H, Dk), std=s, device=device).to(dt)
    k = _normal(gen, (B, T, H, Dk), std=s, device=device).to(dt)
    v = _normal(gen, (B, T, HV, Dv), device=device).to(dt)
    g = _uniform(gen, (B, T, HV, Dk), g_min, 0.0, device=device).to(dt)
    beta = _uniform(gen, (B, T, HV), 0.0, 1.0, device=device).to(dt)
    S0 = (_normal(gen, (B, HV, Dk, Dv), std=w.s0_std, device=device)
          if w.s0_std is not None else None)
    return {"q": q, "k": k, "v": v, "g": g, "beta": beta, "A_log": None,
            "dt_bias": None, "S0": S0}


def decode_state(w: Workload, seed: Optional[int] = None, device="cpu"):
    """Resident fp32 state S [B,HV,Dk,Dv] ~ N(0, s0_std) for a decode workload."""
    gen = torch.Generator(device=device)
    gen.manual_seed((w.seed if seed is None else seed) * 1000003 + 17)
    return _normal(gen, (w.B, w.HV, w.Dk, w.Dv), std=w.s0_std or 0.0, device=device)


def decode_step_inputs(w: Workload, step: int, seed: Optional[int] = None, device="cpu"):
    """Raw inputs of decode step ``step``: q,k [B,H,Dk], v [B,HV,Dv],
    z [B,HV,Dk], beta-logit [B,HV] in w's dtype; A_log [HV] = 0; dt_bias None."""
    gen = torch.Generator(device=device)
    gen.manual_seed((w.seed if seed is None else seed) * 1000003 + 101 + step)
    dt = w.torch_dtype
    B, H, HV, Dk, Dv = w.B, w.H, w.HV, w.Dk, w.Dv
    q = _normal(gen, (B, H, Dk), device=device).to(dt)
    k = _normal(gen, (B, H, Dk), device=device).to(dt)
    v = _normal(gen, (B, HV, Dv), device=device).to(dt)
    z = _normal(gen, (B, HV, Dk), device=device).to(dt)
    beta = _normal(gen, (B, HV), device=device).to(dt)
    A_log = torch.zeros(HV, dtype=torch.float32, device=device)
    return {"q": q, "k": k, "v": v, "g": z, "beta": beta, "A_log": A_log, "dt_bias": None}
